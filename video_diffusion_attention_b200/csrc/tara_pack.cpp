// tara_pack.cpp -- host packer of the per-token metadata of a packed joint sequence.
//
// A shot is packed as an ordered list of segments (text, native Pictures, the output video,
// the selected motion video, audio, other video references).  Video segments are latent frames
// of patches; every patch token of frame f carries the frame's time on the shared 24 fps clock
// ("TARA: Native Temporal Alignment for MiniMax H3 References", "Wiring it": 24 fps on both
// sides; the guide's temporal RoPE origin is aligned to the output clock, so both videos use
// one clock).  Target tokens carry the binding mask weight ("BFS H3 Reference Attention
// Binding (Experimental)", "Inputs you'll set": no mask, one static mask, or one mask per
// prepared shot frame).
#include <cmath>
#include <cstdint>

#include "tara_attn.h"

namespace {

int check_segment(const tara_segment& s) {
  if (s.kind < 0 || s.kind > TARA_SEG_OTHER_VIDEO) return TARA_ERR_SEGMENT;
  if (s.frames < 1 || s.tokens_per_frame < 1) return TARA_ERR_SEGMENT;
  if (s.kind == TARA_SEG_PICTURE && (s.pic < 1 || s.pic > 9)) return TARA_ERR_SEGMENT;
  if (!std::isfinite(s.t0_s) || !std::isfinite(s.frame_dt_s)) return TARA_ERR_SEGMENT;
  const int64_t len = (int64_t)s.frames * s.tokens_per_frame;
  if (s.mask_len < 0) return TARA_ERR_SEGMENT;
  if (s.mask_len != 0) {
    if (s.kind != TARA_SEG_TARGET || s.mask == nullptr) return TARA_ERR_SEGMENT;
    if (s.mask_len != s.tokens_per_frame && s.mask_len != len) return TARA_ERR_SEGMENT;
  }
  return TARA_OK;
}

}  // namespace

extern "C" {

int64_t tara_packed_length(const tara_segment* segs, int32_t n_segs) {
  if (n_segs < 0) return TARA_ERR_SEGMENT;
  if (n_segs > 0 && segs == nullptr) return TARA_ERR_NULL;
  int64_t total = 0;
  for (int32_t i = 0; i < n_segs; ++i) {
    const int rc = check_segment(segs[i]);
    if (rc != TARA_OK) return rc;
    total += (int64_t)segs[i].frames * segs[i].tokens_per_frame;
    if (total > 0x7fffffffLL) return TARA_ERR_TOO_LARGE;
  }
  return total;
}

int tara_pack_token_meta(const tara_segment* segs, int32_t n_segs, uint8_t* seg, float* time_s,
                         uint8_t* pic, float* m, int32_t N) {
  if (!seg || !time_s || !pic || !m) return TARA_ERR_NULL;
  const int64_t total = tara_packed_length(segs, n_segs);
  if (total < 0) return (int)total;
  if (total != (int64_t)N) return TARA_ERR_CAPACITY;
  int64_t k = 0;
  for (int32_t i = 0; i < n_segs; ++i) {
    const tara_segment& s = segs[i];
    const bool target = s.kind == TARA_SEG_TARGET;
    for (int32_t f = 0; f < s.frames; ++f) {
      const float t = (float)(s.t0_s + (double)f * s.frame_dt_s);
      for (int32_t p = 0; p < s.tokens_per_frame; ++p, ++k) {
        seg[k] = (uint8_t)s.kind;
        time_s[k] = t;
        pic[k] = s.kind == TARA_SEG_PICTURE ? (uint8_t)s.pic : 0;
        float w = 1.0f;
        if (target && s.mask_len != 0)
          w = s.mask_len == s.tokens_per_frame ? s.mask[p]
                                               : s.mask[(int64_t)f * s.tokens_per_frame + p];
        m[k] = w;
      }
    }
  }
  return TARA_OK;
}

}  // extern "C"
