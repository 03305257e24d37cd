"""TARA-biased joint self-attention forward for B200 (sm_100a).

The computation (one joint self-attention layer of a reference-to-video diffusion
transformer): plain scaled dot-product attention over the packed joint token sequence, except
that output-video queries attending to the selected motion video's keys lose
min(strength*(max(dt-window,0)/falloff)^2, cap) on the logit ("TARA: Native Temporal
Alignment for MiniMax H3 References", "The temporal rule"), and output-video queries attending
to Picture i gain m*ln(gain_i) ("BFS H3 Reference Attention Binding (Experimental)",
"The exact rule").  Returns O and the per-row log-sum-exp.

All compute runs in libtara_attn.so (C ABI in include/tara_attn.h); this package only
marshals arguments.  Build the library with `python -m video_diffusion_attention_b200.build`.
"""
from ._binding import (  # noqa: F401
    DeviceMeta, HostMeta, TaraError, attn_forward, attn_forward_host, default_params, device_status, load_library,
    make_params, pack_token_meta, packed_length, params_from, prepare_target_mask,
    quantize_qk_int8, selftest_wait, set_kernel_events, SEG_AUDIO, SEG_GUIDE,
    SEG_OTHER_VIDEO, SEG_PICTURE, SEG_TARGET, SEG_TEXT, TARA_BF16, TARA_FP16, TARA_FP32,
)
