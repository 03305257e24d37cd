"""The C ABI from C (no GPU): a small C99 program includes include/tara_attn.h, links
libtara_attn.so and calls the host-only entry points -- defaults, status names, the packer and
the argument checks of the forward -- so the header is valid C and the boundary works without
Python in between."""
import os
import subprocess

import pytest

from video_diffusion_attention_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <math.h>
#include <stdio.h>
#include <string.h>
#include "tara_attn.h"

static int fail(const char* what) { printf("FAIL %s\n", what); return 1; }

int main(void) {
  tara_params p;
  tara_default_params(&p);
  if (p.window != 0.20f || p.falloff != 0.25f || p.strength != 2.0f || p.cap != 6.0f)
    return fail("defaults");
  if (p.n_extra_bindings != 0 || p.qk_int8 != 0 || p.softmax_scale != 0.0f) return fail("defaults2");
  if (strcmp(tara_status_string(TARA_OK), "ok") != 0) return fail("status");

  /* text 3, Picture 2 x 4, target 2 frames x 3 with a static mask, guide 2 x 3 */
  const float mask[3] = {0.25f, 0.5f, 1.0f};
  tara_segment segs[4];
  memset(segs, 0, sizeof(segs));
  segs[0].kind = TARA_SEG_TEXT;    segs[0].frames = 1; segs[0].tokens_per_frame = 3;
  segs[1].kind = TARA_SEG_PICTURE; segs[1].frames = 1; segs[1].tokens_per_frame = 4; segs[1].pic = 2;
  segs[2].kind = TARA_SEG_TARGET;  segs[2].frames = 2; segs[2].tokens_per_frame = 3;
  segs[2].frame_dt_s = 4.0 / 24.0; segs[2].mask = mask; segs[2].mask_len = 3;
  segs[3].kind = TARA_SEG_GUIDE;   segs[3].frames = 2; segs[3].tokens_per_frame = 3;
  segs[3].t0_s = 1.0 / 24.0; segs[3].frame_dt_s = 4.0 / 24.0;
  const int64_t n = tara_packed_length(segs, 4);
  if (n != 19) return fail("length");
  uint8_t seg[19], pic[19];
  float t[19], m[19];
  if (tara_pack_token_meta(segs, 4, seg, t, pic, m, 19) != TARA_OK) return fail("pack");
  if (seg[0] != TARA_SEG_TEXT || seg[3] != TARA_SEG_PICTURE || pic[3] != 2 || pic[0] != 0)
    return fail("roles");
  if (seg[7] != TARA_SEG_TARGET || m[7] != 0.25f || m[11] != 0.5f || m[12] != 1.0f || m[13] != 1.0f)
    return fail("mask");
  if (t[10] != (float)(4.0 / 24.0) || t[13] != (float)(1.0 / 24.0) ||
      t[16] != (float)(1.0 / 24.0 + 4.0 / 24.0))
    return fail("times");
  if (tara_pack_token_meta(segs, 4, seg, t, pic, m, 18) != TARA_ERR_CAPACITY) return fail("capacity");
  segs[1].pic = 10;
  if (tara_packed_length(segs, 4) != TARA_ERR_SEGMENT) return fail("segment");

  /* the forward rejects bad arguments before touching any device */
  if (tara_attn_forward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) != TARA_ERR_NULL)
    return fail("null");
  tara_tensor q = {(void*)0x10000, TARA_BF16, 1, 2, 19, 96};
  tara_token_meta meta;
  memset(&meta, 0, sizeof(meta));
  meta.seg = seg; meta.time_s = t; meta.pic = pic; meta.m = m; meta.N = 19;
  if (tara_attn_forward(&q, &q, &q, &meta, &p, &q, (float*)0x20000, NULL) != TARA_ERR_HEAD_DIM)
    return fail("head dim");
  p.falloff = 0.0f;
  q.D = 128;
  if (tara_attn_forward(&q, &q, &q, &meta, &p, &q, (float*)0x20000, NULL) != TARA_ERR_PARAM)
    return fail("param");
  printf("OK\n");
  return 0;
}
"""


def test_c_program_uses_the_abi(tmp_path):
    lib = libbuild.build()
    src = tmp_path / "caller.c"
    exe = tmp_path / "caller"
    src.write_text(PROGRAM)
    libdir = os.path.dirname(lib)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(exe), "-L", libdir, "-ltara_attn",
                           "-Wl,-rpath," + libdir, "-lm"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "OK", out.stdout + out.stderr
